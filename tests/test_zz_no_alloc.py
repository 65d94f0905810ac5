"""he_rescale_noalloc: the rescale for callers that must not allocate device
memory while they run.  It must give the same residues as he_rescale (the
bit-exact bar of every parity test here), on two calls in a row that share
its fixed scratch array, and must not change the device's free memory: not
on its first call on a freshly created context either (the context's
creation loads its kernels and looks up its array, which CUDA would
otherwise do lazily on first use).

This file is collected last so that a failure here does not stop the rest of
the GPU suite; it also passes when run alone in a fresh process."""
import numpy as np
import pytest
import torch

from oracle import ckks as C
import seeded_inputs as S
from tests.helpers import Setup, lib

pytestmark = pytest.mark.gpu


def _random_ct(P, level, seed):
    c = S.uniform_residues(seed, "ct_residues", P.q[:level], P.N, lead=(2,))
    return C.make_ct(c, level, 2.0 ** 80)


@pytest.mark.parametrize("log_n,L,K,level", [(16, 24, 8, 24), (12, 3, 1, 3), (11, 7, 3, 5)])
def test_noalloc_rescale_matches_he_rescale_twice(log_n, L, K, level):
    he = lib()
    st = Setup(log_n, L, K, 3, seed=900 + log_n)
    P = st.P
    outs = []
    for call in range(2):
        ct = _random_ct(P, level, 1000 * log_n + call)
        x = st.to_gpu(ct)
        y = st.empty_gpu(level)
        # call 0 is the context's first call of any entry point that launches work
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        he.he_rescale_noalloc(st.ctx, x, y)
        he.he_sync(st.ctx)
        assert torch.cuda.mem_get_info()[0] == free_before, call
        ref = st.to_gpu(ct)
        he.he_rescale(st.ctx, ref)  # the existing entry point, in place
        he.he_sync(st.ctx)
        assert y.level == level - 1 and y.scale == ref.scale
        got, want = st.from_gpu(y), st.from_gpu(ref)
        assert np.array_equal(got, want)
        # and the oracle agrees
        assert np.array_equal(got, C.rescale(ct, P)["c"])
        outs.append(got)
    assert not np.array_equal(outs[0], outs[1])


def test_noalloc_rescale_rejects_bad_calls():
    he = lib()
    st = Setup(12, 3, 1, 3, seed=5)
    P = st.P
    x = st.to_gpu(_random_ct(P, 3, 1))
    with pytest.raises(he.HEError) as ei:
        he.he_rescale_noalloc(st.ctx, x, x)  # output overlaps input
    assert ei.value.code == he.HE_EINVAL
    one = st.to_gpu(_random_ct(P, 1, 2))
    y = st.empty_gpu(3)
    with pytest.raises(he.HEError) as ei:
        he.he_rescale_noalloc(st.ctx, one, y)
    assert ei.value.code == he.HE_ELEVEL
