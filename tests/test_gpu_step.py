"""A whole decode step (block install, both views over every layer, consensus,
commit) through the device-resident driver, eager and replayed from CUDA
graphs, against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from lossless_diffusion_speculative_b200 import binding as ob
from lossless_diffusion_speculative_b200 import workloads as wl
from lossless_diffusion_speculative_b200.step import DecodeStep
from gpu_util import assert_attn_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("order,chunk", [("cold", 0), ("interleaved", 0), ("cold", 2), ("cold", (1, 2)),
                                         ("cold", {"diff": (1, 2), "ar": 3})])
@pytest.mark.parametrize("graph", [False, True])
def test_step_matches_oracle(order, chunk, graph):
    # chunk: each view as layer groups (install, then attention, per group),
    # the segmentation the end-to-end benchmark feeds from the host (a group
    # size, or group sizes with the last repeated)
    w = wl.WORKLOADS["qwen3_8b_step"].with_(ctx_lo=1500, ctx_hi=1500, layers=3,
                                            plant="fixed:9")
    st = DecodeStep(w, order=order)
    if graph:
        s = torch.cuda.Stream()
        graphs = st.capture(s, chunk=chunk)
        with torch.cuda.stream(s):
            for _, g in graphs:
                g.replay()
    else:
        st.run_eager(chunk)
    res = st.result()
    assert int(st.status.item()) == 0
    ci = st.consensus_in
    np.testing.assert_array_equal(res.accepted, ci.planted_accept)
    np.testing.assert_array_equal(res.next_token, ci.planted_next)
    np.testing.assert_array_equal(res.ctx_after, w.ctx_lens() + np.minimum(ci.planted_accept + 1, w.K))
    # the last layer's outputs of both views (block of each view installed)
    last = w.layers - 1
    for view in (ob.DIFF, ob.AR):
        li = wl.layer_inputs(w, last, view, poison=False)
        ref = oracle.attention(view, li.q, li.k_cache, li.v_cache, li.ctx_lens)
        assert_attn_close(st.out[view].cpu().numpy(), ref, f"step/{order}/{view}")
