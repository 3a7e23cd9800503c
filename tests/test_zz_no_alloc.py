"""gsq_uniforms_noalloc: the step's Philox uniforms for callers that cannot
call cudaMalloc (their device memory is reserved by another allocator, or
their framework forbids device allocation on its execution path).  Its device
staging is a fixed array inside the library instead of an allocation; this
checks, through the C ABI, that two calls in a row return exactly what the
allocating entry point gsq_debug_uniforms returns (uniforms are bit-exact),
that they equal the oracle's Philox uniforms directly (including counters
whose low word wraps past 2^32), and that counts above the array's capacity
are refused."""
import ctypes as C

import numpy as np
import pytest

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


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_noalloc_uniforms_match_allocating_entry_point(g, mode):
    import torch
    from post_weight_quantization_philox_b200 import synth
    seed = 0x0123_4567_89AB_CDEF
    cfg = synth.small_config(8, 128, 8, mode)
    lay = g.gsq_init(torch.from_numpy(synth.make_weight(cfg)).cuda(),
                     torch.from_numpy(synth.make_calib(cfg)).cuda(), 128, mode,
                     seed=seed)
    L = g.NUM_LOGITS[mode]
    lib = g.lib()
    # two calls in a row; the second is smaller, so stale scratch contents
    # from the first would show up if they leaked into the output
    for t, c0, n in [(3, 1000, g.GSQ_NOALLOC_MAX_COORDS), (9, (1 << 32) - 5, 777)]:
        ref = lay.uniforms(t, c0, n)
        out = np.full((n, L), -1.0, np.float32)
        st = lib.gsq_uniforms_noalloc(mode, seed, t, c0, n, out.ctypes.data, None)
        assert st == g.GSQ_OK, g.error_string(st)
        assert np.array_equal(out.view(np.uint32), ref.view(np.uint32))
    # directly against the oracle's uniforms (the oracle is test
    # infrastructure: plain C from the published Philox definition), across
    # the 2^32 boundary of the counter's low word
    import oracle
    for t, c0, n in [(0, 0, 4096), (12, (1 << 32) - 2048, 4096)]:
        out = np.full((n, L), -1.0, np.float32)
        st = lib.gsq_uniforms_noalloc(mode, seed, t, c0, n, out.ctypes.data, None)
        assert st == g.GSQ_OK, g.error_string(st)
        ref = oracle.uniforms(mode, seed, t, c0, n)
        assert np.array_equal(out.view(np.uint32), ref.view(np.uint32))
    # device output buffer
    dev = torch.zeros((513, L), dtype=torch.float32, device="cuda")
    st = lib.gsq_uniforms_noalloc(mode, seed, 4, 77, 513, dev.data_ptr(), None)
    assert st == g.GSQ_OK
    assert np.array_equal(dev.cpu().numpy().view(np.uint32),
                          lay.uniforms(4, 77, 513).view(np.uint32))
    lay.close()


def test_noalloc_rejects_counts_beyond_capacity(g):
    lib = g.lib()
    out = np.zeros((2, 5), np.float32)
    big = g.GSQ_NOALLOC_MAX_COORDS + 1
    assert lib.gsq_uniforms_noalloc(2, 0, 0, 0, big, out.ctypes.data, None) == g.GSQ_ERR_INVALID_ARG
    assert lib.gsq_uniforms_noalloc(7, 0, 0, 0, 2, out.ctypes.data, None) == g.GSQ_ERR_INVALID_ARG
    assert lib.gsq_uniforms_noalloc(0, 0, 0, 0, 0, out.ctypes.data, None) == g.GSQ_ERR_INVALID_ARG
    assert lib.gsq_uniforms_noalloc(0, 0, 0, 0, 2, None, None) == g.GSQ_ERR_INVALID_ARG
