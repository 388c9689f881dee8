"""Host-side sampler entry points of the C ABI (no GPU needed): the logit-normal
schedule and the guidance schedule against the oracle, and argument checks."""

import numpy as np
import pytest

from oracle import ig4_sampler as S
from tests.gpu_common import lib


@pytest.fixture(scope="module")
def ig4():
    return lib()


@pytest.mark.parametrize("n,mu,std,h,w", [(48, 0.0, 1.5, 1024, 1024), (20, 0.0, 1.75, 512, 512),
                                          (12, 0.5, 1.75, 2048, 352), (1, 0.0, 1.0, 512, 512),
                                          (1000, 0.1, 1.2, 1024, 768), (5, 3.0, 0.3, 256, 256)])
def test_flow_schedule_matches_oracle(ig4, n, mu, std, h, w):
    got = np.array(ig4.ig4_flow_schedule(n, mu, std, h, w))
    ref = S.flow_schedule(n, mu, std, h, w)
    assert got[0] == 1.0 and got[-1] == 0.0
    assert np.max(np.abs(got - ref)) <= 1e-13


@pytest.mark.parametrize("name", sorted(S.PRESETS))
def test_guidance_schedule_presets(ig4, name):
    p = S.PRESETS[name]
    got = ig4.ig4_guidance_schedule(p["num_steps"], p["n_polish"], S.GW_MAIN, S.GW_POLISH)
    assert got == list(S.guidance_schedule(p["num_steps"], p["n_polish"]))


def test_schedule_argument_errors(ig4):
    for args in [(0, 0.0, 1.0, 512, 512), (4, 0.0, 0.0, 512, 512), (4, 0.0, -1.0, 512, 512),
                 (4, float("nan"), 1.0, 512, 512), (4, 0.0, 1.0, 0, 512)]:
        with pytest.raises(ig4.Ig4Error) as e:
            ig4.ig4_flow_schedule(*args)
        assert e.value.status == ig4.IG4_ERR_INVALID_ARG
    with pytest.raises(ig4.Ig4Error) as e:
        ig4.ig4_guidance_schedule(4, 5)
    assert e.value.status == ig4.IG4_ERR_INVALID_ARG
