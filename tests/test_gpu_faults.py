"""Failure handling through the C ABI, without faulting, trapping or hanging
the GPU.

* Allocation failure: the library's pool is told (host side) to fail the
  k-th next allocation, for every k until an init needs fewer; each init
  must return GSQ_ERR_OOM with *out NULL and leave the pool's handed-out
  bytes exactly where they were (nothing leaks on any error path), and a
  clean init must follow.
* Bounded device waits: a context's next forward GEMM is told to wait, with a
  short bound, on a barrier that nothing arrives at, before it issues any
  load or MMA.  The wait runs out; the step must surface GSQ_ERR_TIMEOUT at
  the next sync, the context must then refuse work (sticky GSQ_ERR_STATE),
  and a fresh context on the same device must run a clean step that equals
  an untouched context's.  Needs a B200."""
import ctypes as C

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


def used(g):
    import torch
    b = C.c_uint64()
    assert g.lib().gsq_debug_pool_used(torch.cuda.current_device(), C.byref(b)) == g.GSQ_OK
    return b.value


def every_allocation_fails_cleanly(g, make, limit=200):
    """Fails allocation k of make() for k = 0, 1, ... until make() succeeds;
    returns the number of allocations make() performs."""
    base = used(g)
    try:
        for k in range(limit):
            g.lib().gsq_debug_fail_alloc(k)
            try:
                obj = make()
            except g.GSQError as e:
                assert e.status == g.GSQ_ERR_OOM, (k, e)
                assert used(g) == base, f"allocation {k}: {used(g) - base} bytes leaked"
                continue
            g.lib().gsq_debug_fail_alloc(-1)
            assert k > 0
            obj.close()
            assert used(g) == base
            return k
        raise AssertionError("make() never succeeded")
    finally:
        g.lib().gsq_debug_fail_alloc(-1)


@pytest.mark.parametrize("mode,state16", [(0, False), (2, False), (1, True)])
def test_layer_init_allocation_failures(g, mode, state16):
    import torch
    cfg = synth.small_config(200, 384, 136, mode, number=95)
    W = torch.from_numpy(synth.make_weight(cfg)).cuda()
    X = torch.from_numpy(synth.make_calib(cfg)).cuda()
    n = every_allocation_fails_cleanly(
        g, lambda: g.gsq_init(W, X, 128, mode, seed=1, state_bf16=state16))
    assert n >= 10  # the context's buffers, its staging, the debug words
    # the hook is off again: a normal init and step
    lay = g.gsq_init(W, X, 128, mode, seed=1, state_bf16=state16)
    lay.run(np.array([1.0, 0.5], np.float32), 1e-3)
    assert np.isfinite(lay.last_loss())
    lay.close()


def test_mlp_stage_init_allocation_failures(g):
    import torch
    Xn, Wg, Wu, Wd = synth.make_mlp_stage(128, 256, 384, seed=5)
    R = np.zeros((128, 256), np.float32)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    args = [dev(a) for a in (Xn, R, Wg, Wu, Wd)]
    n = every_allocation_fails_cleanly(g, lambda: g.gsq_mlp_init(*args, grid_mode=0, seed=2))
    assert n >= 10


def test_gptq_workspace_allocation_failure(g):
    import torch
    cfg = synth.small_config(128, 256, 128, 0, number=96)
    W = torch.from_numpy(synth.make_weight(cfg)).cuda()
    X = torch.from_numpy(synth.make_calib(cfg)).cuda()
    base = used(g)
    g.lib().gsq_debug_fail_alloc(0)
    try:
        with pytest.raises(g.GSQError) as e:
            g.gsq_gptq(W, X, 128, 0)
        assert e.value.status == g.GSQ_ERR_OOM
    finally:
        g.lib().gsq_debug_fail_alloc(-1)
    assert used(g) == base
    lev, sc = g.gsq_gptq(W, X, 128, 0)
    assert lev.shape == (128, 256)


def test_bounded_wait_timeout_is_reported_and_sticky(g):
    import torch
    cfg = synth.small_config(256, 512, 256, 0, number=97)
    W = torch.from_numpy(synth.make_weight(cfg)).cuda()
    X = torch.from_numpy(synth.make_calib(cfg)).cuda()
    taus = np.array([1.0, 0.7, 0.5], np.float32)
    ref = g.gsq_init(W, X, 128, 0, seed=4)
    ref.run(taus, 1e-3)
    ref_loss = ref.last_loss()
    ref_logits = ref.get(g.GSQ_DBG_LOGITS)
    ref.close()

    lay = g.gsq_init(W, X, 128, 0, seed=4)
    lay.run(taus[:1], 1e-3)
    assert np.isfinite(lay.last_loss())
    lib = g.lib()
    assert lib.gsq_debug_stall_probe(lay.ctx) == g.GSQ_OK
    # the step itself only enqueues work
    assert lib.gsq_step(lay.ctx, 0.7, 1e-3, 0.9, 0.99) == g.GSQ_OK
    loss = C.c_double()
    assert lib.gsq_last_loss(lay.ctx, C.byref(loss)) == g.GSQ_ERR_TIMEOUT
    # sticky: every later call refuses
    assert lib.gsq_step(lay.ctx, 0.5, 1e-3, 0.9, 0.99) == g.GSQ_ERR_STATE
    assert lib.gsq_last_loss(lay.ctx, C.byref(loss)) == g.GSQ_ERR_STATE
    assert lib.gsq_debug_stall_probe(lay.ctx) == g.GSQ_ERR_STATE
    lay.close()

    # the device is fine: a fresh context follows the untouched one exactly
    again = g.gsq_init(W, X, 128, 0, seed=4)
    again.run(taus, 1e-3)
    assert again.last_loss() == ref_loss
    assert np.array_equal(again.get(g.GSQ_DBG_LOGITS), ref_logits)
    again.close()
