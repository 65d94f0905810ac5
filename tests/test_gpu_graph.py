"""CUDA graph capture of a launch-bound sequence (the tiny configuration,
N = 2^12: NTT round trip, three rotations, one HMult-relin-rescale): the
calls captured on the context's stream and replayed give the eager calls'
residues, and a replay after the input is overwritten in place gives the
oracle's result for the new input.  A call that would grow its scratch
during a capture is refused before any CUDA work."""
import numpy as np
import pytest
import torch

from oracle import ckks as C
import seeded_inputs as S
from tests.helpers import Setup, lib

pytestmark = pytest.mark.gpu

STEPS = (1, 2, -1)


def _sequence(he, ctx, x, d, outs):
    he.he_ntt_inv(ctx, d, 1, 3, 0)
    he.he_ntt_fwd(ctx, d, 1, 3, 0)
    for s_, y in zip(STEPS, outs[:3]):
        he.he_rotate(ctx, x, s_, y)
    he.he_hmult_relin_rescale(ctx, x, x, outs[3])


def test_graph_replay_matches_eager_and_oracle():
    he = lib()
    st = Setup(12, 3, 1, 3, seed=S.master_seed(0))
    P = st.P
    for s_ in STEPS:
        st.upload_rot(s_)
    st.upload_relin()
    z = S.complex_slots(st.seed, P.n_slots, -1, 1)
    ct = st.encrypt(z, 3)
    x = st.to_gpu(ct)
    d = torch.from_numpy(S.uniform_residues(st.seed, "ntt_residues", P.q[:3], P.N).view(np.int64).copy()).cuda()
    d0 = d.clone()

    eager = [st.empty_gpu(3) for _ in range(4)]
    _sequence(he, st.ctx, x, d, eager)  # also sizes the scratch
    he.he_sync(st.ctx)
    assert torch.equal(d, d0)  # NTT round trip

    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    outs = [st.empty_gpu(3) for _ in range(4)]
    g = torch.cuda.CUDAGraph()
    he.he_set_stream(st.ctx, cap)
    with torch.cuda.stream(cap):
        g.capture_begin()
        _sequence(he, st.ctx, x, d, outs)
        g.capture_end()
    he.he_set_stream(st.ctx, torch.cuda.current_stream())
    torch.cuda.current_stream().wait_stream(cap)

    g.replay()
    torch.cuda.synchronize()
    for a, b in zip(outs, eager):
        assert a.level == b.level and a.scale == b.scale
        assert torch.equal(a.data, b.data)
    assert torch.equal(d, d0)

    # a new input written in place: the replay reads it
    z2 = S.complex_slots(st.seed, P.n_slots, -1, 1, 7)
    ct2 = st.encrypt(z2, 3, ct_id=7)
    x.data.copy_(st.to_gpu(ct2).data)
    g.replay()
    torch.cuda.synchronize()
    for s_, y in zip(STEPS, outs[:3]):
        assert np.array_equal(st.from_gpu(y), C.rotate(ct2, s_, st.oracle_rot_key(s_), P)["c"])
    want = C.hmult_relin_rescale(ct2, ct2, st.oracle_relin_key(), P)
    assert np.array_equal(st.from_gpu(outs[3]), want["c"])
    del g


@pytest.mark.filterwarnings("ignore:The CUDA Graph is empty")
def test_capture_refuses_scratch_growth():
    he = lib()
    st = Setup(12, 3, 1, 3, seed=S.master_seed(0))
    st.upload_rot(1)
    x = st.to_gpu(st.encrypt(S.complex_slots(st.seed, st.P.n_slots, -1, 1), 3))
    y = st.empty_gpu(3)
    he.he_sync(st.ctx)
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    he.he_set_stream(st.ctx, cap)
    with torch.cuda.stream(cap):
        g.capture_begin()
        with pytest.raises(he.HEError) as ei:  # no eager run yet: the rotation's scratch would grow
            he.he_rotate(st.ctx, x, 1, y)
        g.capture_end()
    he.he_set_stream(st.ctx, torch.cuda.current_stream())
    assert ei.value.code == he.HE_EINVAL
    assert "capture" in he.he_last_error(st.ctx)
    # outside the capture the same call runs
    he.he_rotate(st.ctx, x, 1, y)
    he.he_sync(st.ctx)
    del g
