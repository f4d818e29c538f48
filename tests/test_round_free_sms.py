"""The round's choice of SMs the draft leaves to the side stream (host logic).

The one-launch draft gives each group of 128 requests (SMs - free) / groups
CTAs, which split the vocabulary's 256-entry tiles; the draft's time follows
the most tiles any CTA streams. The round leaves the most SMs free (up to its
cap) that keep that maximum within 8/7 of the maximum at the library's default
of 2 free SMs."""
import pytest

from speculative_decoding_draft_sample_b200 import spec_round as sr
from speculative_decoding_draft_sample_b200 import workloads as wl


def _brute_tiles(num_sms, B, V, free):
    # every CTA's share, enumerated: CTA c of a group takes tiles c, c + per_m, ...
    m = -(-B // 128)
    n = -(-V // 256)
    free = min(max(free, 0), num_sms - m)
    per_m = max(1, (num_sms - free) // m)
    return max(len(range(c, n, per_m)) for c in range(per_m))


@pytest.mark.parametrize("B,V", [(256, 129280), (64, 151936), (128, 151936), (1024, 151936),
                                 (300, 76760), (4, 1024), (129, 300)])
def test_tiles_per_cta_matches_enumeration(B, V):
    for free in (0, 2, 12, 20, 40, 146, 10000):
        assert sr.draft_tiles_per_cta(148, B, V, free) == _brute_tiles(148, B, V, free), (B, V, free)


def test_choices_at_the_benchmark_shapes():
    # DSpark-5: 505 tiles per group of 128 requests, 73 CTAs per group -> 7 tiles;
    # 20 free SMs -> 64 CTAs -> 8 tiles (8 <= 7 * 8/7)
    assert sr.draft_tiles_per_cta(148, 256, 129280, 2) == 7
    assert sr.beside_free_sms(148, 256, 129280) == 20
    assert sr.draft_tiles_per_cta(148, 256, 129280, 20) == 8
    # one group over V = 151936 (594 tiles): 5 tiles per CTA with 2 or with 29 free
    # (119 CTAs), 6 with 30 free (118 CTAs)
    for B in (64, 128):
        assert sr.beside_free_sms(148, B, 151936) == 29
        assert sr.draft_tiles_per_cta(148, B, 151936, 29) == 5
        assert sr.draft_tiles_per_cta(148, B, 151936, 30) == 6
    # Stress: 8 groups, 18 CTAs each -> 33 tiles; 12 free -> 17 CTAs -> 35 <= 37;
    # 13 free -> 16 CTAs -> 38 > 37
    assert sr.beside_free_sms(148, 1024, 151936) == 12
    assert sr.draft_tiles_per_cta(148, 1024, 151936, 13) == 38


@pytest.mark.parametrize("w", list(wl.ALL.values()), ids=lambda w: w.name)
def test_choice_is_within_the_slack_and_the_cap(w):
    f = sr.beside_free_sms(148, w.B, w.V)
    assert sr.DEFAULT_FREE_SMS <= f <= sr.MAX_FREE_SMS
    t0 = sr.draft_tiles_per_cta(148, w.B, w.V, sr.DEFAULT_FREE_SMS)
    assert sr.draft_tiles_per_cta(148, w.B, w.V, f) <= t0 * sr.FREE_SMS_SLACK + 1e-9
    # no larger count within the cap keeps the bound
    for g in range(f + 1, sr.MAX_FREE_SMS + 1):
        assert sr.draft_tiles_per_cta(148, w.B, w.V, g) > t0 * sr.FREE_SMS_SLACK + 1e-9
