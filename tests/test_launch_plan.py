"""The sampler's launch planning on the host (no device): which scheme a batch
gets, the cluster sizes and parts of both kernels, and the grid of the pass
over marked rows, through ``vsl_sample_plan_for``."""
import pytest

import vocab_sharded_logits_b200 as vsl

PREFERRED_PART, MAX_PART = 20480, 32768


def _expected(R, V, sms, maxc):
    c = 1
    while c < 16 and -(-V // c) > PREFERRED_PART:
        c *= 2
    while c > maxc:
        c //= 2
    part = -(-(-(-V // c)) // 4) * 4
    sc = max([x for x in (1, 2, 4, 8) if R * x <= 2 * sms] or [1])
    side = R <= sms
    return {
        "launches": 3 if side else 2, "side_by_side": int(side),
        "stream_cluster": sc, "stream_part": -(-(-(-V // sc)) // 4) * 4, "stream_grid": R * sc,
        "cluster": c, "part": part, "others_grid": R * c if side else 0,
        "deferred_grid": max(1, min(R, 2 * sms // c)) * c,
    }


@pytest.mark.parametrize("R", [1, 8, 64, 74, 148, 149, 512, 9600])
@pytest.mark.parametrize("S,V_s", [(4, 37984), (8, 31040), (8, 32768), (8, 18992), (2, 512)])
@pytest.mark.parametrize("sms,maxc", [(148, 16), (148, 8), (132, 8)])
def test_plan_matches_the_rules(R, S, V_s, sms, maxc):
    V = S * V_s
    got = vsl.sample_plan(R, S, V_s, sms, maxc)
    assert got == _expected(R, V, sms, maxc)
    # what the rules are for
    assert got["cluster"] * got["part"] >= V and got["part"] % 4 == 0 and got["part"] <= MAX_PART
    assert got["stream_cluster"] * got["stream_part"] >= V
    assert got["deferred_grid"] <= max(2 * sms, got["cluster"])
    if got["side_by_side"]:
        assert got["stream_cluster"] >= 2 and got["stream_grid"] <= 2 * sms
    else:
        assert got["stream_cluster"] == 1  # one CTA per row: the streaming kernel also takes top-k-off rows


def test_the_configurations_on_a_148_sm_part():
    decode = vsl.sample_plan(64, 4, 37984, 148, 16)
    assert decode["launches"] == 3 and decode["stream_cluster"] == 4 and decode["cluster"] == 8
    assert decode["part"] == 18992 and decode["deferred_grid"] == 296
    spec = vsl.sample_plan(512, 4, 37984, 148, 16)
    assert spec["launches"] == 2 and spec["stream_grid"] == 512 and spec["deferred_grid"] == 296
    wide = vsl.sample_plan(64, 8, 31040, 148, 16)
    assert wide["cluster"] == 16 and wide["part"] == 15520 and wide["deferred_grid"] == 18 * 16
    assert vsl.sample_plan(64, 8, 31040, 148, 8)["part"] == 31040


@pytest.mark.parametrize("args,status", [
    ((0, 4, 1024, 148, 8), "VSL_ERR_INVALID_ARG"),
    ((4, 0, 1024, 148, 8), "VSL_ERR_INVALID_ARG"),
    ((4, 4, 1024, 0, 8), "VSL_ERR_INVALID_ARG"),
    ((4, 4, 1024, 148, 0), "VSL_ERR_INVALID_ARG"),
    ((4, 4, 1022, 148, 8), "VSL_ERR_ALIGNMENT"),
    ((4, 17, 1024, 148, 8), "VSL_ERR_UNSUPPORTED"),
    ((4, 16, 65536, 148, 16), "VSL_ERR_UNSUPPORTED"),   # 2^20 logits: more than 16 parts of 32,768
    ((4, 16, 32768, 148, 8), "VSL_ERR_UNSUPPORTED"),    # 2^19 logits on clusters of at most 8
])
def test_plan_rejects_what_vsl_sample_rejects(args, status):
    with pytest.raises(vsl.VslError) as e:
        vsl.sample_plan(*args)
    assert status in str(e.value)
