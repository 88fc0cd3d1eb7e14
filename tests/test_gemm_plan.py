"""owq_gemm_plan, the prefill product's launch shape, on the host (no GPU needed).

The plan is a model, so these tests pin what holds for any sensible choice -- token tile
widths, every split non-empty with at least 4 steps, no tail when the last wave of whole tiles
is (nearly) full, a tail where it is short -- plus the choices on the LLaMA-13B layer pair that
bench.py times."""
import itertools

import pytest

from tests.test_abi import owq  # noqa: F401  (module fixture: builds and loads the library)

SMS = 148   # B200


def _plan(owq, N, K, M, sms=SMS):
    st, p = owq.owq_gemm_plan(N, K, M, sms)
    assert st == 0, (N, K, M, sms)
    return p


def test_errors(owq):
    assert owq.owq_gemm_plan(0, 128, 1, SMS)[0] == 2          # N < 1
    assert owq.owq_gemm_plan(128, 100, 1, SMS)[0] == 2        # K not a multiple of 128
    assert owq.owq_gemm_plan(128, 65536 + 128, 1, SMS)[0] == 2
    assert owq.owq_gemm_plan(128, 128, 0, SMS)[0] == 2        # M < 1
    assert owq.owq_gemm_plan(128, 128, 65537, SMS)[0] == 2
    assert owq.owq_gemm_plan(128, 128, 1, 0)[0] == 12         # sms < 1
    assert owq.LIB.owq_gemm_plan(128, 128, 1, SMS, None) == 1  # OWQ_ERR_NULL


def test_tile_width(owq):
    for M, bn in ((1, 64), (64, 64), (65, 128), (256, 128), (257, 256), (65536, 256)):
        assert _plan(owq, 4096, 4096, M)["tile_tokens"] == bn


@pytest.mark.parametrize("N,K", [(128, 128), (4096, 4096), (5120, 13824), (13824, 5120), (2816, 4096),
                                 (5100, 4096), (131072, 128), (40, 65536)])
def test_invariants(owq, N, K):
    nK = K // 128
    for M, sms in itertools.product((1, 17, 64, 100, 256, 300, 1000, 2048, 4096, 65536), (1, 16, 132, 148)):
        p = _plan(owq, N, K, M, sms)
        bn = p["tile_tokens"]
        tiles = -(-N // 128) * -(-M // bn)
        assert p["splits"] == 1 or p["tail_tiles"] == 0    # never both
        if tiles >= sms:
            assert p["splits"] == 1
        for sp in (p["splits"], p["tail_splits"]):
            assert 1 <= sp <= max(1, nK // 4)
            if sp > 1:                                      # the splits formed, each at least 4 steps
                ks = -(-nK // sp)
                assert -(-nK // ks) == sp and ks >= 4
        if p["tail_tiles"]:
            assert p["tail_splits"] > 1 and tiles > sms
            assert 1 <= p["tail_tiles"] < -(-M // bn)
            assert tiles % sms != 0                         # whole waves leave nothing idle
        else:
            assert p["tail_splits"] == 1


def test_few_tiles_split_every_tile(owq):
    p = _plan(owq, 5120, 13824, 64)        # 40 tiles on 148 SMs
    assert p["splits"] == 3 and p["tail_tiles"] == 0
    p = _plan(owq, 128, 128, 1)            # one step of K: nothing to split
    assert p["splits"] == 1


def test_tail_where_the_last_wave_is_short(owq):
    # LLaMA-13B down 5120 x 13824 at 2048 tokens: 40 x 8 = 320 tiles = 2 waves + 24 tiles
    p = _plan(owq, 5120, 13824, 2048)
    assert p["tail_tiles"] == 1 and p["tail_splits"] >= 2
    # LLaMA-13B up 13824 x 5120: 864 tiles = 5 waves + 124 (the last wave 84% full): unsplit
    p = _plan(owq, 13824, 5120, 2048)
    assert p["tail_tiles"] == 0 and p["splits"] == 1
    # exact waves: 148 x 2 tiles
    p = _plan(owq, 148 * 128, 4096, 512)
    assert p["tail_tiles"] == 0
