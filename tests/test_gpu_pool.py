"""The library's device memory pool (gsq_pool.cu): contexts built in memory
that an earlier context freed, or after the reserve went back to the driver,
behave exactly like the first one.  Needs a B200."""
import numpy as np
import pytest

from post_weight_quantization_philox_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from post_weight_quantization_philox_b200 import build
    build.build()
    from post_weight_quantization_philox_b200 import gsq
    return gsq


def trajectory(g, W, X, mode, taus):
    import torch
    lay = g.gsq_init(torch.from_numpy(W).cuda(), torch.from_numpy(X).cuda(), 128, mode, seed=7)
    lay.run(taus, 1e-3)
    out = [lay.get(w) for w in (g.GSQ_DBG_LOGITS, g.GSQ_DBG_MOM, g.GSQ_DBG_SCALES)]
    out.append(lay.last_loss())
    return lay, out


@pytest.mark.parametrize("mode", [0, 2])
def test_reused_and_released_memory(g, mode):
    cfg = synth.small_config(256, 512, 192, mode, number=95, outlier_cols=4, outlier_scale=10.0)
    W, X = synth.make_weight(cfg), synth.make_calib(cfg)
    taus = synth.tau_schedule(1.0, 0.05, 8)
    a, ra = trajectory(g, W, X, mode, taus)
    # a second context while the first is alive, then one in the first's memory
    b, rb = trajectory(g, W, X, mode, taus)
    a.close()
    c, rc = trajectory(g, W, X, mode, taus)
    b.close()
    c.close()
    g.gsq_release_cached_memory()
    d, rd = trajectory(g, W, X, mode, taus)
    d.close()
    # with no reserve kept, every context maps fresh memory
    g.gsq_set_cached_memory_limit(0)
    try:
        e, re_ = trajectory(g, W, X, mode, taus)
        e.close()
        f, rf = trajectory(g, W, X, mode, taus)
        f.close()
    finally:
        g.gsq_set_cached_memory_limit(2 ** 64 - 1)
    for other in (rb, rc, rd, re_, rf):
        for x, y in zip(ra, other):
            assert np.array_equal(np.asarray(x), np.asarray(y))
