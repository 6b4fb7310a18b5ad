"""The allocation-free timestep entry point (h3dit_time_embed_static) gives the
same result as the context-based one (h3dit_time_embed).

Some callers cannot allocate device memory at all (a plugin that may only touch
the buffers its host application hands it, or a serving process that forbids
allocation after start-up), so they cannot lend a context its workspace; this
entry point keeps its scratch in a fixed array inside the library instead. The
test calls it twice in a row through the C ABI, each time against the
workspace-based entry point on the same inputs, and checks that sizes past the
array are refused before anything runs. It passes on its own in a fresh
process as well as after the other tests.
"""
import ctypes as C

import pytest

from image_generation_b200 import synth
from oracle import dit_block as O
from tests.helpers import assert_close, time_tensors, to_np

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.mark.parametrize("dims", [synth.SMALL, synth.FULL_96], ids=["hidden768", "hidden5376"])
def test_static_time_embed_matches_context_entry_point(dims):
    from image_generation_b200 import h3dit as H

    tw_np = synth.time_weights(dims, 21)
    tw = time_tensors(tw_np)
    bw = {k: torch.zeros(16, device="cuda", dtype=torch.bfloat16) for k in
          ("w_qkv", "w_o", "w_ff1", "w_ff2", "w_ada")}
    bw["b_ada"] = torch.zeros(16, device="cuda")
    cfg = H.make_config(dims.hidden, dims.heads, dims.head_dim, dims.ffn, 1, 16)
    ctx = H.Context(cfg, tw, [bw])
    stream = torch.cuda.current_stream().cuda_stream
    D = dims.hidden
    for t in (0.25, 0.8):  # two calls in a row on the shared scratch array
        want = torch.empty(D, device="cuda")
        got = torch.full((D,), float("nan"), device="cuda")
        ctx.time_embed(t, want)
        st = H.lib.h3dit_time_embed_static(tw["w_t1"].data_ptr(), tw["b_t1"].data_ptr(),
                                           tw["w_t2"].data_ptr(), tw["b_t2"].data_ptr(), D, t,
                                           cfg.t_scale, got.data_ptr(), stream)
        assert st == H.H3DIT_OK
        torch.cuda.synchronize()
        assert ctx.sync_status() == 0
        assert_close(to_np(got), to_np(want), f"static vs context time embed, t={t}",
                     cos_min=0.999999, rel_max=1e-4)
        ocfg = O.config_for(D, dims.heads, dims.head_dim, dims.ffn)
        assert_close(to_np(got), O.timestep_condition(t, tw_np, ocfg), "static time embed vs oracle",
                     cos_min=0.999999, rel_max=1e-4)
    ctx.close()


def test_static_time_embed_refuses_sizes_past_its_scratch():
    from image_generation_b200 import h3dit as H

    big = H.H3DIT_STATIC_TIME_MAX_HIDDEN
    buf = torch.zeros(64, device="cuda")
    p = buf.data_ptr()
    stream = torch.cuda.current_stream().cuda_stream
    assert H.lib.h3dit_time_embed_static(p, p, p, p, big + 4, 0.5, 1000.0, p, stream) \
        == H.H3DIT_ERR_UNSUPPORTED
    assert H.lib.h3dit_time_embed_static(p, p, p, p, 6, 0.5, 1000.0, p, stream) \
        == H.H3DIT_ERR_INVALID_ARG
    assert H.lib.h3dit_time_embed_static(None, p, p, p, 64, 0.5, 1000.0, p, stream) \
        == H.H3DIT_ERR_INVALID_ARG
    torch.cuda.synchronize()
